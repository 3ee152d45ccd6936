import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: oracle-heavy CPU work (full-size parity)")


def read_golden(name):
    """Parse a `key = value` fixture; '#' starts a comment."""
    out = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line or "=" not in line:
                continue
            k, v = line.split("=", 1)
            out[k.strip()] = v.strip()
    return out


def floats(s):
    return [float(t) for t in s.replace(";", " ").split()]


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


def cuda_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def qlib():
    """The CUDA library through its Python binding; GPU tests only."""
    if not cuda_available():
        pytest.skip("no CUDA device")
    import bit_nf4_quantized_22_b200 as q
    q.load()
    return q
