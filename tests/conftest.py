import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size checks (minutes)")


def dense_mask_eventwise(events, b, N):
    """Visibility written straight from the replay rule, one event at a time:
    start from the causal mask and, for every event of sequence b, hide its
    range from every query at or after its time. Independent of the oracle's
    kill-time formulation."""
    m = np.tril(np.ones((N, N), dtype=bool))
    for (s, tau, a, e) in np.asarray(events).reshape(-1, 4):
        if s == b:
            m[tau:, a:e] = False
    return m


def pytest_terminal_summary(terminalreporter):
    """Parity report of the GPU comparisons: per check family the largest flat
    max |got - want| next to the largest excess beyond the stored value's
    rounding (what the assertions bound). Also written as JSON lines to
    $KVS_PARITY_REPORT when that is set."""
    gu = sys.modules.get("gpu_util")
    if gu is None or not gu.REPORT:
        return
    fam = {}
    for what, flat, exc, tol in gu.REPORT:
        # one row per check family and tolerance (bf16 and fp32 runs of a check apart)
        key = (what.split(" b")[0].split(" call")[0], tol)
        f0, e0, n0 = fam.get(key, (0.0, -1e30, 0))
        fam[key] = (max(f0, flat), max(e0, exc), n0 + 1)
    tr = terminalreporter
    tr.write_sep("-", "parity: flat max-abs | excess beyond rounding | tolerance (checks)")
    for key in sorted(fam):
        f, e, n = fam[key]
        tr.write_line(f"{key[0][:48]:48s} {f:10.3g} {e:10.3g} {key[1]:8.2g} ({n})")
    path = os.environ.get("KVS_PARITY_REPORT")
    if path:
        import json
        with open(path, "w") as fh:
            for what, flat, exc, tol in gu.REPORT:
                fh.write(json.dumps({"check": what, "flat_max_abs": flat, "excess": exc, "tol": tol}) + "\n")


@pytest.fixture
def rng():
    return np.random.default_rng(1234)
