"""Shared pytest configuration: the ``gpu`` marker and common helpers."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an NVIDIA B200 (sm_100a) GPU")


def golden_path(name: str) -> str:
    return os.path.join(ROOT, "tests", "golden", name)


def read_golden_numbers(name: str):
    vals = []
    with open(golden_path(name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                vals.extend(line.split())
    return vals


@pytest.fixture(scope="session")
def gpu_lib():
    """The CUDA library, built in-tree; fails loudly when it is missing."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_fully_quantized_b200 as F
    F.load()
    return F
