import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def build_lib():
    """Builds libspx.so in-tree (without importing the package, which needs it)."""
    import importlib.util
    path = os.path.join(ROOT, "long_context_decode_indexpool_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_spx_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session")
def golden_constants():
    path = os.path.join(ROOT, "tests", "golden", "page_constants.txt")
    out = {}
    with open(path, encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs = line.split("|", 1)[0]
            k, v = lhs.split("=")
            out[k.strip()] = int(v.strip())
    return out
