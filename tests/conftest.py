import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")
    config.addinivalue_line("markers", "slow: CPU test that takes more than a few seconds")


@pytest.fixture(scope="session")
def toy():
    import gen
    return gen.workload_inputs("toy")


def _numpy_oracle():
    """The numpy oracle under the names the C++ oracle's wrapper uses."""
    from types import SimpleNamespace
    from oracle import e4m3, moe
    ns = SimpleNamespace(**{k: getattr(moe, k) for k in dir(moe) if not k.startswith("_")})
    ns.e4m3_table = lambda: e4m3.DECODE
    ns.e4m3_decode = e4m3.decode
    ns.e4m3_encode = e4m3.encode
    ns.name = "numpy"
    return ns


def _cpp_oracle():
    from oracle import cpp
    cpp.name = "cpp"
    return cpp


@pytest.fixture(scope="session", params=["numpy", "cpp"])
def O(request):
    """Each oracle pin runs on both oracle implementations: the numpy one and
    the plain-loop C++ one."""
    return _numpy_oracle() if request.param == "numpy" else _cpp_oracle()
