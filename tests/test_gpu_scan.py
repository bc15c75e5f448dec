"""GPU parity of the chunked SSD scan (and of the full prefill layer) against
the fp64 oracle on identical seeded inputs, called through the C ABI.

Sizes span several chunks and a ragged last chunk; the full-size workloads
are checked element by element (configs 0-2) or on a 4096-token prefix plus
size-independent properties (the 262144-token one).  Both tensor-core
kernels are covered: dense batches whose groups hold an even number of
heads run head pairs (e.g. 2, 4, 6, 8 and 16 heads per group below, the
8B and long-context workloads), the others one head per item (1, 3 and 5
heads per group, the 3B workload); each in its dense and long-chain forms,
with long-memory heads (|A| down to 0.01) and with strong decay (|A| up to
50, dt up to 2.1), where the decay factors of masked-out columns overflow."""
import math

import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_output, assert_state, cuda, f64, norm_max_abs
from ssd_selective_scan_b200 import layer, synth

pytestmark = pytest.mark.gpu


def _oracle_scan(inp, s, L=None):
    L = s.L if L is None else L
    x, B, C = synth.split_channels(inp["u"][:, :L], s)
    return oracle.selective_scan(
        f64(x).reshape(s.b, L, s.H, s.P), f64(B).reshape(s.b, L, s.G, s.N),
        f64(C).reshape(s.b, L, s.G, s.N), f64(inp["dt_raw"][:, :L]), f64(inp["A"]),
        f64(inp["dt_bias"]), f64(inp["D"]),
        None if inp["init_state"] is None else f64(inp["init_state"]))


def _gpu_scan(inp, s, u=None, L=None, init_state="inp", final_state=True):
    L = s.L if L is None else L
    # the ABI takes one token stride and batch stride L * row_stride
    ud = cuda(inp["u"][:, :L]) if u is None else u.contiguous()
    x, B, C = layer.split_channels(ud, s.H, s.P, s.G, s.N)
    init = cuda(inp["init_state"]) if isinstance(init_state, str) else init_state
    dt = cuda(inp["dt_raw"][:, :L].contiguous())
    y, fs = layer.chunk_scan_fwd(x, B, C, dt, cuda(inp["A"]), cuda(inp["dt_bias"]),
                                 cuda(inp["D"]), init, Q=s.Q, final_state=final_state)
    return y, fs


def _check(y, fs, y_ref, fs_ref, s, what):
    torch.cuda.synchronize()
    e = assert_output(y, y_ref, s.dtype, f"{what} y")
    es = assert_state(fs, fs_ref, s.dtype, f"{what} final state")
    return e, es


CASES = {
    "tiny_fp32": (synth.CONFIGS[0], {}),
    "f32_ragged_n128": (synth.CONFIGS[0].with_(b=2, L=200, H=4, N=128, G=2), dict(init_state=True)),
    "bf16_ragged_q128": (synth.CONFIGS[1].with_(b=2, L=300, H=8, G=2), dict(init_state=True)),
    "bf16_q64_g_eq_h": (synth.CONFIGS[1].with_(b=1, L=200, H=4, G=4, Q=64), {}),
    # the tensor-core path (bf16, P 64, N 128, Q 128) with one head per group
    # and with two: every head runs its own recurrence on its group's B and C
    "bf16_tc_g_eq_h": (synth.CONFIGS[1].with_(b=2, L=300, H=8, G=8), dict(init_state=True)),
    "bf16_tc_two_heads_per_group": (synth.CONFIGS[1].with_(b=2, L=300, H=8, G=4), dict(dt_bias=True)),
    "bf16_g1": (synth.CONFIGS[1].with_(b=1, L=256, H=6, G=1), dict(dt_bias=True)),
    "bf16_long_memory": (synth.CONFIGS[1].with_(b=1, L=640, H=4, G=2),
                         dict(a_range=(0.01, 2.0), init_state=True)),
    "bf16_short_L": (synth.CONFIGS[1].with_(b=3, L=5, H=4, G=2), dict(init_state=True)),
    "bf16_n16": (synth.CONFIGS[1].with_(b=1, L=130, H=4, N=16, G=1), {}),
    # more (sequence, head) chains than the persistent grid has CTAs: chains
    # are cut between CTAs and finished from a handed-over state
    "bf16_many_chains_handoff": (synth.CONFIGS[1].with_(b=3, L=300, H=128, G=8), dict(init_state=True)),
    "bf16_many_chains_long_memory": (synth.CONFIGS[1].with_(b=5, L=520, H=64, G=8),
                                     dict(a_range=(0.01, 2.0))),
    # strong decay (|A| 12 to 50, dt 0.7 to 2.1: the state keeps between
    # 2^-12 and 2^-153 of itself per token), so the decay factors of
    # masked-out columns overflow and those of early columns underflow; head
    # pairs and one head per item
    "bf16_tc_strong_decay_pairs": (synth.CONFIGS[1].with_(b=2, L=300, H=8, G=4),
                                   dict(a_range=(8.0, 64.0), dt_range=(0.0, 2.0), init_state=True)),
    "bf16_tc_strong_decay_one_head": (synth.CONFIGS[1].with_(b=2, L=300, H=6, G=2),
                                      dict(a_range=(8.0, 64.0), dt_range=(0.0, 2.0), init_state=True)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_scan_matches_oracle(name):
    s, kw = CASES[name]
    inp = synth.scan_inputs(s, 31000 + len(name), **kw)
    y_ref, fs_ref = _oracle_scan(inp, s)
    y, fs = _gpu_scan(inp, s)
    _check(y, fs, y_ref, fs_ref, s, name)


@pytest.mark.parametrize("cfg", [0, 1, 2])
def test_scan_full_size_matches_oracle(cfg):
    s = synth.CONFIGS[cfg]
    inp = synth.scan_inputs(s, synth.config_seed(cfg))
    y_ref, fs_ref = _oracle_scan(inp, s)
    y, fs = _gpu_scan(inp, s)
    _check(y, fs, y_ref, fs_ref, s, s.name)


def test_long_context_prefix_causality_and_handoff():
    """262144 tokens: the oracle checks a 4096-token prefix (y and state from a
    separate 4096-token call); the full call must reproduce that prefix's y
    bit for bit (causality, same chunking: no range of the full call starts
    inside its first 4096 tokens), two sampled heads of the full call match
    the oracle over all 262144 tokens (the full call cuts every chain into
    ranges that rebuild their starting states), and a hand-off at token
    131072 through init_state must reproduce the full call's second half."""
    s = synth.CONFIGS[3]
    inp = synth.scan_inputs(s, synth.config_seed(3))
    Lp = 4096
    y_ref, fs_ref = _oracle_scan(inp, s, L=Lp)
    ud = cuda(inp["u"])
    yp, fsp = _gpu_scan(inp, s, u=ud[:, :Lp], L=Lp)
    _check(yp, fsp, y_ref, fs_ref, s.with_(L=Lp), "prefix")
    y, fs = _gpu_scan(inp, s, u=ud)
    torch.cuda.synchronize()
    assert torch.equal(y[:, :Lp], yp), "full call's prefix differs from the prefix call"
    # heads 5 and 42 (groups 0 and 5) over the whole sequence, one by one
    heads, hpg = [5, 42], s.H // s.G
    x, B, C = synth.split_channels(inp["u"], s)
    x = x.reshape(s.b, s.L, s.H, s.P)[:, :, heads]
    B = B.reshape(s.b, s.L, s.G, s.N)[:, :, [h // hpg for h in heads]]
    C = C.reshape(s.b, s.L, s.G, s.N)[:, :, [h // hpg for h in heads]]
    ys_ref, fss_ref = oracle.selective_scan(
        f64(x), f64(B), f64(C), f64(inp["dt_raw"][:, :, heads]), f64(inp["A"][heads]),
        f64(inp["dt_bias"][heads]), f64(inp["D"][heads]), None)
    del x, B, C
    _check(y[:, :, heads], fs[:, heads], ys_ref, fss_ref, s, "sampled heads, full length")
    half = s.L // 2
    _, f_half = _gpu_scan(inp, s, u=ud[:, :half], L=half)
    inp2 = dict(inp, dt_raw=inp["dt_raw"][:, half:])
    y2, fs2 = _gpu_scan(inp2, s.with_(L=s.L - half), u=ud[:, half:], init_state=f_half)
    torch.cuda.synchronize()
    assert norm_max_abs(y2, y[:, half:]) <= 1e-2
    assert norm_max_abs(fs2, fs) <= 1e-3
    assert torch.isfinite(y).all()


LONG = {
    # fewer chains than SMs: each chain is cut into equal ranges of >= 32
    # chunks, and each range after the first rebuilds its starting state
    # from the 32 chunks before it (2 chains of 157 chunks -> 4 ranges each)
    "rebuilt_start": (synth.CONFIGS[1].with_(b=1, L=20000, H=2, G=1), dict(init_state=True)),
    # 2 chains of 64 chunks -> 2 ranges each: the second starts at chunk 32,
    # so its walk back reaches the chain's start and adds the decayed
    # initial state
    "walk_reaches_chain_start": (synth.CONFIGS[1].with_(b=1, L=8100, H=2, G=2),
                                 dict(init_state=True, dt_bias=True)),
    # long-memory heads (|A| down to 0.01): over 32 chunks their decay stays
    # above 2^-64, so those ranges wait for the state published before them;
    # the other heads rebuild theirs
    "long_memory_falls_back": (synth.CONFIGS[1].with_(b=2, L=30000, H=4, G=2),
                               dict(a_range=(0.01, 2.0), init_state=True)),
    # 32 chains of 256 chunks (32 heads in 4 groups): 4 aligned ranges per
    # chain, 128 CTAs, with an initial state and dt_bias
    "aligned_ranges_32_heads": (synth.CONFIGS[1].with_(b=1, L=32768, H=32, G=4),
                                dict(init_state=True, dt_bias=True)),
    # head pairs (2 heads per group): 2 pair chains of 64 chunks -> 2 ranges
    # each; the second range's walk reaches the chain's start and adds both
    # heads' decayed initial states
    "pairs_walk_reaches_chain_start": (synth.CONFIGS[1].with_(b=1, L=8100, H=4, G=2),
                                       dict(init_state=True, dt_bias=True)),
    # one head per item (3 heads per group) with long-memory heads: 6 chains
    # of 157 chunks, 4 ranges each, some rebuilt and some waiting for the
    # published state
    "odd_groups_long_memory": (synth.CONFIGS[1].with_(b=1, L=20000, H=6, G=2),
                               dict(a_range=(0.01, 2.0), init_state=True)),
    # head pairs with strong decay: every rebuilding walk stops after its
    # first chunk, whose decay already falls below 2^-64 for both heads
    "pairs_strong_decay_cut": (synth.CONFIGS[1].with_(b=1, L=8100, H=4, G=2),
                               dict(a_range=(8.0, 64.0), dt_range=(0.0, 2.0), init_state=True)),
}


@pytest.mark.parametrize("name", sorted(LONG))
def test_long_chains_match_oracle(name):
    s, kw = LONG[name]
    inp = synth.scan_inputs(s, 61000 + len(name), **kw)
    y_ref, fs_ref = _oracle_scan(inp, s)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ud = cuda(inp["u"])
    x, B, C = layer.split_channels(ud, s.H, s.P, s.G, s.N)
    y, fs = layer.chunk_scan_fwd(x, B, C, cuda(inp["dt_raw"]), cuda(inp["A"]), cuda(inp["dt_bias"]),
                                 cuda(inp["D"]), cuda(inp["init_state"]), Q=s.Q, status=status)
    _check(y, fs, y_ref, fs_ref, s, name)
    assert int(status.item()) == 0, "a bounded wait gave up"


def test_split_prefill_and_decode_extend_prefill():
    """prefill(0..t) then prefill(t..L) from its state, and prefill(L-1) then a
    decode step, agree with one prefill(L) and with the oracle."""
    s = synth.CONFIGS[1].with_(b=2, L=385, H=8, G=2)
    inp = synth.scan_inputs(s, 555, init_state=True)
    y_ref, fs_ref = _oracle_scan(inp, s)
    ud = cuda(inp["u"])
    t = 200
    ya, fa = _gpu_scan(inp, s.with_(L=t), u=ud[:, :t], L=t)
    inp_b = dict(inp, dt_raw=inp["dt_raw"][:, t:])
    yb, fb = _gpu_scan(inp_b, s.with_(L=s.L - t), u=ud[:, t:], init_state=fa)
    _check(torch.cat([ya, yb], 1), fb, y_ref, fs_ref, s, "split prefill")
    L1 = s.L - 1
    _, f1 = _gpu_scan(inp, s.with_(L=L1), u=ud[:, :L1], L=L1)
    xd, Bd, Cd = layer.split_channels(ud[:, L1], s.H, s.P, s.G, s.N)
    yd = layer.state_update(f1, xd, Bd, Cd, cuda(inp["dt_raw"][:, L1].contiguous()),
                            cuda(inp["A"]), cuda(inp["dt_bias"]), cuda(inp["D"]))
    torch.cuda.synchronize()
    assert norm_max_abs(yd, y_ref[:, L1]) <= 2e-2
    assert norm_max_abs(f1, fs_ref) <= 2e-2


def test_empty_sequence_copies_state():
    s = synth.CONFIGS[1].with_(b=2, L=0, H=8, G=2)
    init = torch.randn(2, 8, 64, 128, device="cuda")
    x = torch.zeros(2, 0, s.conv_dim, dtype=torch.bfloat16, device="cuda")
    xv, Bv, Cv = layer.split_channels(x, s.H, s.P, s.G, s.N)
    dt = torch.zeros(2, 0, 8, dtype=torch.bfloat16, device="cuda")
    A = -torch.ones(8, device="cuda")
    y, fs = layer.chunk_scan_fwd(xv, Bv, Cv, dt, A, init_state=init)
    torch.cuda.synchronize()
    assert y.numel() == 0 and torch.equal(fs, init)


def test_layer_prefill_matches_oracle():
    """conv1d+SiLU then the scan, against the oracle run from the raw xBC
    (so the bf16 rounding of the conv output is inside the bound too)."""
    s = synth.CONFIGS[1].with_(b=2, L=520)
    inp = synth.layer_inputs(s, 777, conv_bias=True, conv_state=True, init_state=True)
    y_ref, fs_ref, cs_ref = oracle.layer_prefill(
        f64(inp["xBC"]), f64(inp["w"]), f64(inp["bias"]), f64(inp["conv_state"]),
        f64(inp["dt_raw"]), f64(inp["A"]), f64(inp["dt_bias"]), f64(inp["D"]),
        f64(inp["init_state"]), s.H, s.P, s.G, s.N)
    cs = cuda(inp["conv_state"])
    y, fs = layer.layer_prefill(cuda(inp["xBC"]), cuda(inp["w"]), cuda(inp["dt_raw"]),
                                cuda(inp["A"]), s.H, s.P, s.G, s.N, bias=cuda(inp["bias"]),
                                conv_state=cs, dt_bias=cuda(inp["dt_bias"]), D=cuda(inp["D"]),
                                init_state=cuda(inp["init_state"]), Q=s.Q)
    _check(y, fs, y_ref, fs_ref, s, "layer prefill")
    assert np.array_equal(f64(cs), cs_ref)


def test_scan_is_deterministic():
    s = synth.CONFIGS[1].with_(b=2, L=512, H=16)
    inp = synth.scan_inputs(s, 99)
    y1, f1 = _gpu_scan(inp, s)
    y2, f2 = _gpu_scan(inp, s)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(f1, f2)
