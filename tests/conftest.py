import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")


_CACHE = {}


@pytest.fixture(scope="session")
def inputs_cache():
    """Session cache of seeded inputs: key (config, experts) -> dict of arrays."""
    import workloads

    def get(cfg, experts=True):
        key = (cfg, experts)
        if key not in _CACHE:
            if (cfg, True) in _CACHE:
                return _CACHE[(cfg, True)]
            _CACHE[key] = workloads.make_inputs(cfg, experts=experts)
        return _CACHE[key]

    return get
