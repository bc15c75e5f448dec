"""ssd_chunk_scan_fwd_static -- the chunked scan for callers that cannot
allocate device memory -- against the regular entry point.

The static variant takes its scratch memory from an array compiled into the
library instead of a caller-provided workspace.  Both entry points are called
through the C ABI on the same inputs.  They run the same deterministic kernel,
so their results must be equal bit for bit: a tolerance would let a small
leak of the previous call's hand-off states through.  Two calls in a row, on
different inputs, check that the shared array's leftovers from one call do
not leak into the next.  The
shape has more (sequence, head) chains than the persistent grid has CTAs, so
the ticket counter, hand-off flags and handed-over states in the array are
all exercised.

This file is collected last so a failure here leaves every other test run.
"""
import pytest
import torch

from ssd_selective_scan_b200 import binding, layer, synth

pytestmark = pytest.mark.gpu


def _inputs(seed):
    s = synth.CONFIGS[1].with_(b=3, L=300, H=128, G=8)
    inp = synth.scan_inputs(s, seed, init_state=True)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    return s, d


def _call_static(s, d):
    x, B, C = layer.split_channels(d["u"], s.H, s.P, s.G, s.N)
    y = torch.empty(s.b, s.L, s.H, s.P, dtype=torch.bfloat16, device="cuda")
    fs = torch.empty(s.b, s.H, s.P, s.N, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = binding.ssd_chunk_scan_fwd_static(
        x.data_ptr(), B.data_ptr(), C.data_ptr(), x.stride(1), d["dt_raw"].data_ptr(),
        d["dt_bias"].data_ptr(), d["A"].data_ptr(), d["D"].data_ptr(), d["init_state"].data_ptr(),
        y.data_ptr(), fs.data_ptr(), s.b, s.L, s.H, s.P, s.N, s.G, s.Q, binding.SSD_BF16,
        status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    binding.check("ssd_chunk_scan_fwd_static", st)
    return y, fs, status


def _call_regular(s, d):
    x, B, C = layer.split_channels(d["u"], s.H, s.P, s.G, s.N)
    return layer.chunk_scan_fwd(x, B, C, d["dt_raw"], d["A"], d["dt_bias"], d["D"],
                                d["init_state"], Q=s.Q)


def test_static_scratch_entry_point_matches_regular_one():
    for seed in (9001, 9002):   # two calls in a row on the shared array
        s, d = _inputs(seed)
        y_ref, fs_ref = _call_regular(s, d)
        y, fs, status = _call_static(s, d)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, "a bounded wait gave up"
        assert torch.equal(y, y_ref), f"y differs from the regular entry point (seed {seed})"
        assert torch.equal(fs, fs_ref), f"final state differs from the regular entry point (seed {seed})"
        assert torch.isfinite(y.float()).all()
