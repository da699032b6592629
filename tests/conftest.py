import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _ensure_built():
    """Build the generator, the oracle and the CUDA library if they are missing or stale."""
    import importlib.util
    import seeded_inputs
    import oracle
    seeded_inputs.build()
    oracle.build()
    spec = importlib.util.spec_from_file_location(
        "na_build", os.path.join(ROOT, "neighborhood_attention_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


_ensure_built()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on CPU")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.load()
