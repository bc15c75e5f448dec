"""Write the oracle regression fixtures in this folder.

Calls only ``oracle`` (and fixed literal inputs), so every stored value comes
from the fp64 oracle, whose arithmetic is pinned by tests/oracle_checks.py.
The fixtures then guard the oracle against silent drift: a later change to its
arithmetic must regenerate them, and its commit must say why.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def tiny_layer_case():
    """One small layer call: conv1d(k=4)+SiLU over x|B|C, then the scan.
    Recurrence: "Hybrid Architectures for Language Models" summary page,
    section 2 Background; conv over x, B and C with a k-column cache: the same
    page, appendix C (Mamba cache size)."""
    rng = np.random.default_rng(20260099)
    b, L, H, P, N, G, k = 1, 9, 2, 2, 3, 1, 4
    cd = H * P + 2 * G * N
    inp = {
        "xBC": np.round(rng.standard_normal((b, L, cd)), 3),
        "w": np.round(rng.standard_normal((cd, k)) * 0.5, 3),
        "bias": np.round(rng.standard_normal(cd) * 0.3, 3),
        "conv_state": np.round(rng.standard_normal((b, cd, k)), 3),
        "dt_raw": np.round(rng.uniform(-4, 1, (b, L, H)), 3),
        "dt_bias": np.round(rng.standard_normal(H) * 0.5, 3),
        "A": np.round(-np.exp(rng.uniform(0, np.log(16), H)), 3),
        "D": np.round(rng.standard_normal(H), 3),
        "init_state": np.round(rng.standard_normal((b, H, P, N)) * 0.3, 3),
    }
    y, fs, cs = oracle.layer_prefill(inp["xBC"], inp["w"], inp["bias"], inp["conv_state"],
                                     inp["dt_raw"], inp["A"], inp["dt_bias"], inp["D"],
                                     inp["init_state"], H, P, G, N, nthreads=1)
    return {
        "citation": tiny_layer_case.__doc__.strip(),
        "shape": dict(b=b, L=L, H=H, P=P, N=N, G=G, k=k),
        "inputs": {k_: v.tolist() for k_, v in inp.items()},
        "expected": {"y": y.tolist(), "final_state": fs.tolist(), "conv_state_out": cs.tolist()},
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_tiny_layer.json"), "w") as f:
        json.dump(tiny_layer_case(), f, indent=1)
    print("wrote oracle_tiny_layer.json")
