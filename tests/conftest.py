import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a B200)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle_mod():
    mutant = os.environ.get("QMM_ORACLE_MUTANT_SRC")
    if mutant:
        # tests/test_oracle_mutations.py: the pins run against a copy of the oracle's C source
        # with one planted mistake, built beside that copy (a separate module instance)
        import importlib.util
        spec = importlib.util.spec_from_file_location("oracle_mutant", os.path.join(ROOT, "oracle", "__init__.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod._SRC = mutant
        mod._LIB_PATH = os.path.splitext(mutant)[0] + ".so"
        mod._lib = None
        mod.build(force=True)
        return mod
    import oracle
    oracle.build()
    return oracle
