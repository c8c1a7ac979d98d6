import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload parity (minutes)")


def ensure_built():
    """Build libsage.so if a source is newer (loads build.py by path, so the
    package, which loads the library, is not imported first)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_sage_build", os.path.join(ROOT, "action_diffusion_transformers_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="session")
def adt():
    """The CUDA library binding; it raises ImportError when libsage.so is missing."""
    ensure_built()
    import action_diffusion_transformers_b200 as m
    return m
