import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: multi-GB layer shapes")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def moe():
    """The CUDA library's binding, for GPU tests (fails when there is no device)."""
    import torch
    import top_routing_grouped_03_b200 as m
    m.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def golden(name: str) -> dict:
    """Parse a ``key = value  # comment`` fixture from tests/golden/."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name), encoding="utf-8") as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line or "=" not in line:
                continue
            k, v = line.split("=", 1)
            out[k.strip()] = v.strip()
    return out


def size_bytes(text: str) -> float:
    num, unit = text.split()
    return float(num) * {"B": 1, "KiB": 2 ** 10, "MiB": 2 ** 20, "GiB": 2 ** 30}[unit]
