import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: longer CPU test")


@pytest.fixture(scope="session")
def oracle():
    import oracle as _oracle
    _oracle.build()
    return _oracle


@pytest.fixture(autouse=True)
def _checks_build_sites(request):
    """Under the checks build (DFW_LIBRARY=checks), every GPU test also fails
    if any range check of the kernels fired while it ran."""
    yield
    if os.environ.get("DFW_LIBRARY", "") != "checks" or request.node.get_closest_marker("gpu") is None:
        return
    import ctypes

    import lossless_entropy_coded_canonical_b200 as dfw
    enabled, site = ctypes.c_uint32(0), ctypes.c_uint32(0)
    assert dfw.lib().dfw_checks_report(ctypes.byref(enabled), ctypes.byref(site)) == dfw.OK
    assert enabled.value == 1, "DFW_LIBRARY=checks but the library has no checks"
    assert site.value == 0, f"a range check failed at site {site.value}"
