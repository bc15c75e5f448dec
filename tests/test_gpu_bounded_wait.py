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

from parity_util import TOL_BF16_NMA, norm_max_abs
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
    y2, _ = layer.chunk_scan_fwd(x, B, C, d["dt_raw"], d["A"], d["dt_bias"], d["D"], None, Q=s.Q)
    assert norm_max_abs(y, y2) <= TOL_BF16_NMA
    assert torch.isfinite(y.float()).all()
