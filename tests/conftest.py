import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: large host-side work (full-size workloads)")


@pytest.fixture(scope="session")
def oracle():
    import oracle as o
    o.lib()
    return o


_PROBLEMS = {}


@pytest.fixture(scope="session")
def problem_cache():
    """Seeded workloads are costly to draw at full size; share them across tests."""
    from synth import make_problem

    def get(name, **kw):
        key = (name, tuple(sorted(kw.items())))
        if key not in _PROBLEMS:
            _PROBLEMS[key] = make_problem(name, **kw)
        return _PROBLEMS[key]
    return get


@pytest.fixture(scope="session")
def qgmm():
    """The binding over the in-tree CUDA library (built here if missing or stale)."""
    from quantized_moe_grouped_persistent_b200 import build
    build.build()
    import quantized_moe_grouped_persistent_b200 as q
    q.lib()
    return q
