"""Failure detection on the GPU without a fault: a bounded wait runs out.

Every device wait of the tensor-core scan gives up after a time limit,
records SSD_ERR_TIMEOUT in the call's status word and lets its kernel run to
the end.  ssd_selftest_bounded_wait makes that wait run out on purpose (a
barrier nothing arrives on, 5 ms limit).  The test checks the reported
status, that the second wait after the give-up did not wait again (the
self-test reports SSD_ERR_CUDA otherwise), and that the context is still
usable: a scan launched right after gives the oracle's result.
"""
import pytest
import torch

import oracle
from parity_util import assert_output, assert_state, f64
from ssd_selective_scan_b200 import binding, layer, synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = binding.ssd_selftest_bounded_wait(status.data_ptr(), 5_000_000,
                                           torch.cuda.current_stream().cuda_stream)
    binding.check("ssd_selftest_bounded_wait", st)
    torch.cuda.synchronize()
    assert int(status.item()) == binding.SSD_ERR_TIMEOUT

    # the same context runs a normal scan afterwards, with a clean status
    s = synth.CONFIGS[1].with_(b=1, L=256, H=8, G=2)
    inp = synth.scan_inputs(s, 77)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    x, B, C = layer.split_channels(d["u"], s.H, s.P, s.G, s.N)
    status.zero_()
    y, fs = layer.chunk_scan_fwd(x, B, C, d["dt_raw"], d["A"], d["dt_bias"], d["D"], None, Q=s.Q,
                                 status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    xo, Bo, Co = synth.split_channels(inp["u"], s)
    y_ref, fs_ref = oracle.selective_scan(
        f64(xo).reshape(s.b, s.L, s.H, s.P), f64(Bo).reshape(s.b, s.L, s.G, s.N),
        f64(Co).reshape(s.b, s.L, s.G, s.N), f64(inp["dt_raw"]), f64(inp["A"]), f64(inp["dt_bias"]),
        f64(inp["D"]), None)
    assert_output(y, y_ref, s.dtype, "scan after the self-test: y")
    assert_state(fs, fs_ref, s.dtype, "scan after the self-test: final state")
