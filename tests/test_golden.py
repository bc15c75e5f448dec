"""Oracle regression fixtures (tests/golden/, written by make_golden.py from
the oracle alone) still reproduce: guards the pinned oracle against drift."""
import json
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_tiny_layer_fixture_reproduces():
    with open(os.path.join(GOLDEN, "oracle_tiny_layer.json")) as f:
        fx = json.load(f)
    s = fx["shape"]
    i = {k: np.asarray(v, dtype=np.float64) for k, v in fx["inputs"].items()}
    y, fs, cs = oracle.layer_prefill(i["xBC"], i["w"], i["bias"], i["conv_state"], i["dt_raw"],
                                     i["A"], i["dt_bias"], i["D"], i["init_state"],
                                     s["H"], s["P"], s["G"], s["N"], nthreads=1)
    e = fx["expected"]
    np.testing.assert_allclose(y, e["y"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(fs, e["final_state"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(cs, e["conv_state_out"], rtol=0, atol=0)
