import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_cases(name):
    """Parse a golden file of 'case', then tagged lines of numbers."""
    cases, cur = [], None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tag, _, rest = line.partition(" ")
            if tag == "case":
                cur = {"name": rest}
                cases.append(cur)
            else:
                cur[tag] = np.array([float(v) for v in rest.split()], dtype=np.float64)
    return cases


@pytest.fixture(scope="session")
def c0_layer():
    """Workload c0 (T=64, d=256, h=128) quantised by the oracle's Eq. (6)."""
    import oracle
    from moe_ffn_layer_fp32_b200 import synth
    w = synth.WORKLOADS["c0"]
    lw = synth.workload_layer(w)
    q = oracle.quantize_layer(lw)
    x = synth.workload_x(w)
    return w, lw, q, x


@pytest.fixture(scope="session")
def c0_oracle(c0_layer):
    import oracle
    w, lw, q, x = c0_layer
    y, dumps = oracle.moe_layer(q, x, dumps=True, partials=True)
    return y, dumps
