import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_sessionstart(session):
    # Build the oracle (gcc) and the CUDA library (nvcc cross-compiles without
    # a GPU) if they are missing or older than their sources.
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_nvfp4_build", os.path.join(ROOT, "nvfp4_block_scaled_21_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import oracle
    oracle.build()


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="session")
def facts(golden_dir):
    """Format facts the pages state (tests/golden/format_facts.json, each with its citation)."""
    import json
    with open(os.path.join(golden_dir, "format_facts.json")) as f:
        return json.load(f)


def has_gpu() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False
