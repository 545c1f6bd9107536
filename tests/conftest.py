import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100) GPU")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle.get()


@pytest.fixture(autouse=True)
def _debug_build_checks(request):
    """Under W4_LIBRARY=debug (the index-checking library), every GPU test
    must leave the device error word clear: a failed device-side index check
    records W4_ERR_BOUNDS there."""
    yield
    if os.environ.get("W4_LIBRARY") != "debug" or request.node.get_closest_marker("gpu") is None:
        return
    from w4_quant_matmul_b200 import _lib
    assert _lib.LIB_PATH.endswith("libw4_debug.so")
    rc = _lib.load().w4_check_device_error()
    assert rc == _lib.W4_OK, _lib.status_string(rc)

