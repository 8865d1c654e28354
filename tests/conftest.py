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


@pytest.fixture
def rng():
    return np.random.default_rng(1234)
