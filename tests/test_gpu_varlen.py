"""Ragged prefill (ssd_chunk_scan_fwd_varlen) on the GPU against the oracle.

Sequences of unequal lengths are packed along the token dimension, each
scanned from its own initial state ("Hybrid Architectures for Language
Models", section 2: every sequence is its own recurrence; the serving
reading is a prefill batch of unequal prompts).  The oracle runs each
sequence alone in fp64 on the exact values the GPU consumed.

Covered: the tensor-core path (bf16, P = 64, N = 128, Q = 128) and the
general path (fp32); empty sequences inside and at the end of the batch;
lengths 1, 127/128/129 around a chunk; strong decay; the benchmark's prompt-length
mix; many short sequences (many chains,
tails of 1 token); one long sequence next to short ones, so that scheduling
ranges start and end inside one chain; equal lengths, which must give the
dense call's result bit for bit where both calls take the one-head kernel
(an odd number of heads per group; with an even number the dense call runs
head pairs, whose y is summed in another order, and the two agree within
the bf16 bound); a prompt prefilled as two calls with the
state handed over; and an invalid cu_seqlens, which must write nothing and
report SSD_ERR_INVALID_ARG.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import TOL_BF16_NMA, assert_output, f64, norm_max_abs
from ssd_selective_scan_b200 import binding, layer, synth

pytestmark = pytest.mark.gpu


def _ragged(shape, lens, seed, init=True, dt_bias=True, **decay):
    """Packed inputs of a ragged batch: x [T, H, P], B, C [T, G, N] (views of
    one [T, conv_dim] tensor), dt_raw [T, H], cu_seqlens, per-sequence init.
    dt_bias ~ N(0, 0.5) exercises the bias; dt_bias=False is the workloads'
    recipe (bias 0), which keeps the fp32 cumulative decays in the range the
    1e-4 bound is set for.  `decay` passes a_range / dt_range on."""
    T = int(sum(lens))
    s = shape.with_(b=1, L=max(T, 1))
    inp = synth.scan_inputs(s, seed, dt_bias=dt_bias, **decay)
    u = inp["u"][0, :T].cuda()
    x = u[:, : s.H * s.P].view(T, s.H, s.P)
    B = u[:, s.H * s.P: s.H * s.P + s.G * s.N].view(T, s.G, s.N)
    C = u[:, s.H * s.P + s.G * s.N:].view(T, s.G, s.N)
    dt = inp["dt_raw"][0, :T].contiguous().cuda()
    g = torch.Generator().manual_seed(seed + 1)
    h0 = (torch.randn(len(lens), s.H, s.P, s.N, generator=g) * 0.3).cuda() if init else None
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    return s, dict(x=x, B=B, C=C, dt_raw=dt, A=inp["A"].cuda(), dt_bias=inp["dt_bias"].cuda(),
                   D=inp["D"].cuda(), init_state=h0, cu=cu)


def _run(s, d, **kw):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y, fs = layer.chunk_scan_fwd_varlen(d["x"], d["B"], d["C"], d["dt_raw"], d["A"], d["cu"], d["dt_bias"], d["D"],
                                        d["init_state"], Q=s.Q, status=status, **kw)
    torch.cuda.synchronize()
    return y, fs, int(status.item())


def _oracle(d):
    return oracle.selective_scan_varlen(f64(d["x"]), f64(d["B"]), f64(d["C"]), f64(d["dt_raw"]), f64(d["A"]),
                                        d["cu"].cpu().numpy(), f64(d["dt_bias"]), f64(d["D"]),
                                        None if d["init_state"] is None else f64(d["init_state"]))


def _check(s, d, y, fs, status, dtype):
    assert status == 0
    y_ref, fs_ref = _oracle(d)
    cu = d["cu"].cpu().numpy()
    for i in range(len(cu) - 1):
        a, b = int(cu[i]), int(cu[i + 1])
        if b > a:
            assert_output(y[a:b], y_ref[a:b], dtype, f"y of sequence {i} (length {b - a})")
        # final states: normalised max-abs, as in the dense parity tests
        tol = 1e-4 if dtype == "f32" else TOL_BF16_NMA
        es = norm_max_abs(fs[i], fs_ref[i])
        assert es <= tol, f"final state of sequence {i}: {es:.3e} > {tol}"


BF16 = synth.CONFIGS[1].with_(H=8, G=2)          # tensor-core path: P 64, N 128, Q 128
F32 = synth.CONFIGS[0].with_(H=4, G=2, N=16)     # general path: fp32, Q 64


def test_varlen_tensor_core_path():
    lens = [300, 1, 128, 0, 129, 513, 127, 0]
    s, d = _ragged(BF16, lens, 501)
    y, fs, st = _run(s, d)
    _check(s, d, y, fs, st, "bf16")


def test_varlen_general_path_f32():
    lens = [100, 0, 1, 64, 65, 200, 0]
    s, d = _ragged(F32, lens, 502, dt_bias=False)
    y, fs, st = _run(s, d)
    _check(s, d, y, fs, st, "f32")


def test_varlen_many_short_sequences():
    rng = np.random.default_rng(503)
    lens = list(rng.integers(0, 8, size=300))
    s, d = _ragged(BF16, lens, 503)
    y, fs, st = _run(s, d)
    _check(s, d, y, fs, st, "bf16")


def test_varlen_strong_decay():
    # |A| 12 to 50 and dt 0.7 to 2.1 (no bias): each token keeps between
    # 2^-12 and 2^-153 of the state, so masked-out decay factors overflow
    # and early columns underflow, in full and partial chunks
    lens = [300, 1, 129, 0, 257]
    s, d = _ragged(BF16, lens, 505, dt_bias=False, a_range=(8.0, 64.0), dt_range=(0.0, 2.0))
    y, fs, st = _run(s, d)
    _check(s, d, y, fs, st, "bf16")


def test_varlen_prompt_length_mix():
    # the benchmark's recipe of prompt lengths (log-uniform 64-4096 tokens)
    lens = synth.ragged_lengths(6000, 77)
    assert len(lens) > 2
    s, d = _ragged(BF16, lens, 506)
    y, fs, st = _run(s, d)
    _check(s, d, y, fs, st, "bf16")


def test_varlen_ranges_inside_one_chain():
    # 2 heads x (157 + 1 + 1) chunks over 9 CTAs (fewer chains than SMs, so
    # the long chains are split): ranges start and end inside one chain and
    # rebuild their starting states from the chunks before them
    lens = [20000, 5, 7]
    s, d = _ragged(BF16.with_(H=2, G=1), lens, 504)
    y, fs, st = _run(s, d)
    _check(s, d, y, fs, st, "bf16")


@pytest.mark.parametrize("hpg", [3, 4], ids=["one_head_kernel", "head_pairs"])
def test_varlen_equal_lengths_match_the_dense_call(hpg):
    b, L = 3, 300
    s, d = _ragged(BF16.with_(H=2 * hpg, G=2), [L] * b, 505)
    y, fs, st = _run(s, d)
    assert st == 0
    yd, fsd = layer.chunk_scan_fwd(d["x"].view(b, L, s.H, s.P), d["B"].view(b, L, s.G, s.N),
                                   d["C"].view(b, L, s.G, s.N), d["dt_raw"].view(b, L, s.H), d["A"],
                                   d["dt_bias"], d["D"], d["init_state"], Q=s.Q)
    torch.cuda.synchronize()
    if hpg % 2:   # the same kernel on both calls
        assert torch.equal(y.view(b, L, s.H, s.P), yd)
        assert torch.equal(fs, fsd)
    else:         # the dense call runs head pairs
        assert norm_max_abs(y.view(b, L, s.H, s.P), yd) <= TOL_BF16_NMA
        assert norm_max_abs(fs, fsd) <= TOL_BF16_NMA


def test_varlen_chunked_prefill_hands_the_state_over():
    L, t = 700, 333
    s, d = _ragged(BF16, [L], 506)
    y, fs, _ = _run(s, d)
    first = dict(d, x=d["x"][:t], B=d["B"][:t], C=d["C"][:t], dt_raw=d["dt_raw"][:t].contiguous(),
                 cu=torch.tensor([0, t], dtype=torch.int32, device="cuda"))
    ya, fa, _ = _run(s, first)
    second = dict(d, x=d["x"][t:], B=d["B"][t:], C=d["C"][t:], dt_raw=d["dt_raw"][t:].contiguous(),
                  cu=torch.tensor([0, L - t], dtype=torch.int32, device="cuda"), init_state=fa)
    yb, fb, _ = _run(s, second)
    assert norm_max_abs(torch.cat([ya, yb]), y) <= TOL_BF16_NMA
    assert norm_max_abs(fb, fs) <= TOL_BF16_NMA


@pytest.mark.parametrize("bad", [[0, 50, 40, 100], [1, 50, 100], [0, 50, 99]], ids=["decreasing", "start", "end"])
def test_varlen_invalid_cu_seqlens_writes_nothing(bad):
    s, d = _ragged(BF16, [50, 50], 507)
    d["cu"] = torch.tensor(bad, dtype=torch.int32, device="cuda")
    nseq = len(bad) - 1
    if nseq != 2:
        d["init_state"] = None
    y = torch.full((100, s.H, s.P), 7.0, dtype=torch.bfloat16, device="cuda")
    fs = torch.full((nseq, s.H, s.P, s.N), 7.0, dtype=torch.float32, device="cuda")
    _, _, st = _run(s, d, y=y, final_state=fs)
    assert st == binding.SSD_ERR_INVALID_ARG
    assert bool((y == 7.0).all()) and bool((fs == 7.0).all())
