import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session")
def orc():
    from oracle import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _checked_build_status(request):
    """Under the bounds-checked debug build (NVFP4_LIB=.../libnvfp4_checked.so) every GPU test must
    leave the binding's own status words at 0: no kernel access outside its buffer was skipped
    (and no data-dependent error went unnoticed in a call made without a status argument)."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import bit_kv_cache_24_b200 as nv
    if nv._lib is None or not nv.checked_build():
        return
    code = nv.checked_status()
    assert code == 0, f"checked build: device status {code} ({nv.lib().nvfp4_status_string(code).decode()})"
