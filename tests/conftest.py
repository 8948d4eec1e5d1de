import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


def pytest_collection_modifyitems(config, items):
    # Files named test_zz_* run last so that a run that stops at the first
    # failure has already executed everything else.
    items.sort(key=lambda it: 1 if os.path.basename(str(it.fspath)).startswith("test_zz_") else 0)


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _debug_bounds_sweep(request):
    """With GDN2_DEBUG_BOUNDS=1 every library call goes through the debug build
    (libgdn2_debug.so, device-side range checks); after each GPU test no check
    may have failed.  `GDN2_DEBUG_BOUNDS=1 pytest -m gpu` sweeps the whole suite."""
    yield
    if os.environ.get("GDN2_DEBUG_BOUNDS") != "1" or request.node.get_closest_marker("gpu") is None:
        return
    import gated_delta_rule_92_b200 as g
    assert os.path.basename(g.lib()._name) == "libgdn2_debug.so"
    site = g.debug_bounds_site()
    assert site is None, f"a device-side range check failed: buffer {site[0]}, line {site[1]}"
