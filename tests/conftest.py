import os
import sys

import pytest

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if REPO not in sys.path:
    sys.path.insert(0, REPO)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def built():
    """Builds libmedusa_b200.so and the generator library in-tree (no-op when fresh)."""
    return load_build_module().build_all()


def load_build_module():
    """The build script, loaded by path (the package itself refuses to import
    until the library it builds exists)."""
    import importlib.util
    path = os.path.join(REPO, "speculative_decoding_heads_b200", "_build.py")
    spec = importlib.util.spec_from_file_location("medusa_b200_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod
